"""Sequence-sharded (context-parallel) attention: a ring of K/V chunks.

"【词汇专栏】FlashAttention：大模型训练的加速器" (section 3.2, item 2) splits a
long sequence across devices, each working on its own part, and joins the
parts' attention results.  Adding those results, as the page puts it, is not
attention; the exact join is the log-sum-exp merge of partial results
(fa_lse_merge in include/fa.h), and that is what is done here.

Layout ("zigzag").  With R ranks the sequence of N rows is cut into 2R equal
chunks of C = N / (2R) rows; rank r holds chunks r and 2R-1-r, stored as one
tensor [2, B, H, C, D] (a "shard", chunk r first).  Under causal masking each
rank then owns the same amount of work: one early and one late chunk.

Forward on rank r.  For s = 0 .. R-1 the rank holds the K/V shard of rank
src = (r - s) mod R.  Each of its query chunks a meets each key chunk b of
that shard: b < a is a full (unmasked) square attention, b == a the causal
diagonal, b > a is skipped (non-causal attention takes every pair).  Every
pair is one fa_fwd_merge call on (C x C) chunks, which folds the pair's
(O, LSE) into the query chunk's running fp32 result in its epilogue.  While step s computes, the shard for step
s+1 is already travelling: each rank sends what it holds to rank r+1 and
receives from rank r-1 (NCCL send/recv over NVLink on GPUs, gloo on CPU).

Backward on rank r.  The same pairs, each against the query chunk's FULL
output and LSE (so every pair's dQ, dK, dV are exact terms of the
whole-sequence gradient): the row statistics of each query chunk are formed
once (fa_bwd_stats), and every pair is one fa_bwd_accumulate call that adds
its dQ into the chunk's local fp32 sum and its dK, dV into the fp32 sums of
the K/V shard it holds.  Those sums travel with the shard around the ring and,
after R hops, reach their owner complete.  The next step's K/V transfer
overlaps the current step's kernels; the incoming dK/dV sums are waited for
before the step's pairs add into them.

The per-pair arithmetic, the merge and the accumulation run in the sm_100a
kernels of the C ABI (KernelOps); this module only plans the pairs and moves
chunks.  ``ops`` can be replaced (the tests drive the same schedule with
float64 reference arithmetic on CPU); there is no fallback when it is not.
"""
from __future__ import annotations

import functools
import math
from typing import Sequence

import torch
import torch.distributed as dist


# ------------------------------------------------------------------ layout
def zigzag_chunk_ids(rank: int, world: int) -> tuple[int, int]:
    """The two sequence chunks (of 2 * world) that `rank` holds, early one first."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank, 2 * world - 1 - rank


def chunk_len(N: int, world: int) -> int:
    if N % (2 * world) != 0:
        raise ValueError(f"sequence length {N} must be a multiple of 2 * world = {2 * world}")
    return N // (2 * world)


def shard_sequence(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """[B, H, N, ...] -> this rank's zigzag shard [2, B, H, C, ...] (contiguous)."""
    C = chunk_len(x.shape[2], world)
    a, b = zigzag_chunk_ids(rank, world)
    return torch.stack([x[:, :, a * C:(a + 1) * C], x[:, :, b * C:(b + 1) * C]]).contiguous()


def unshard_sequence(shards: Sequence[torch.Tensor]) -> torch.Tensor:
    """Inverse of shard_sequence over all ranks' shards, in rank order."""
    world = len(shards)
    pieces = [None] * (2 * world)
    for r, s in enumerate(shards):
        a, b = zigzag_chunk_ids(r, world)
        pieces[a], pieces[b] = s[0], s[1]
    return torch.cat(pieces, dim=2)


def pair_plan(rank: int, src: int, world: int, causal: bool) -> list[tuple[int, int, bool]]:
    """(query slot, key slot, causal flag) of every chunk pair that rank `rank`
    computes while it holds the K/V shard of rank `src`; slots index the
    shards' first dimension."""
    qa = zigzag_chunk_ids(rank, world)
    kb = zigzag_chunk_ids(src, world)
    plan = []
    for qs in (0, 1):
        for ks in (0, 1):
            a, b = qa[qs], kb[ks]
            if not causal:
                plan.append((qs, ks, False))
            elif b < a:
                plan.append((qs, ks, False))
            elif b == a:
                plan.append((qs, ks, True))
    return plan


def ring_plans(rank: int, world: int, causal: bool) -> list[tuple[int, list[tuple[int, int, bool]]]]:
    """[(src, pairs)] for steps s = 0 .. world-1 of rank `rank`."""
    out = []
    for s in range(world):
        src = (rank - s) % world
        out.append((src, pair_plan(rank, src, world, causal)))
    return out


def pair_flops(C: int, D: int, B: int, Hq: int, causal_flag: bool, backward: bool) -> float:
    """Flops of one chunk pair under the usual convention: 4 C^2 D per head
    forward, 10 C^2 D backward, half on the causal diagonal."""
    f = (10.0 if backward else 4.0) * C * C * D * B * Hq
    return f / 2 if causal_flag else f


# ------------------------------------------------------------------ arithmetic
class KernelOps:
    """Per-pair arithmetic through the C ABI's sm_100a kernels."""

    acc_dtype = torch.float32

    def __init__(self):
        from . import attention as A  # loads libfa_sm100.so; raises when it is missing
        self.A = A
        self._ws = None

    def empty_acc(self, shape, like: torch.Tensor) -> torch.Tensor:
        return torch.empty(shape, dtype=self.acc_dtype, device=like.device)

    def fwd(self, q, k, v, causal_flag: bool, scale: float):
        return self.A.fwd(q, k, v, causal=causal_flag, scale=scale)

    def bwd(self, q, k, v, o, do, lse, causal_flag: bool, scale: float):
        B, Hq, N, D = q.shape
        need = self.A.workspace_bytes(B, Hq, k.shape[1], N, D, causal_flag, scale)
        if self._ws is None or self._ws.numel() < need or self._ws.device != q.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        return self.A.bwd(q, k, v, o, do, lse, causal=causal_flag, scale=scale, workspace=self._ws)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first: bool, out=None):
        self.A.lse_merge(o_acc, lse_acc, o_part, lse_part, first=first, out=out)

    def fwd_merge(self, q, k, v, causal_flag: bool, scale: float, o_acc, lse_acc, first: bool, out=None):
        self.A.fwd_merge(q, k, v, o_acc, lse_acc, causal=causal_flag, scale=scale, first=first, out=out)

    def bwd_prepare(self, o, do, lse, scale: float):
        return self.A.bwd_stats(o, do, lse, scale=scale)

    def bwd_accumulate(self, q, k, v, do, prep, causal_flag: bool, scale: float, dq_acc, dk_acc, dv_acc,
                       first_dq: bool, first_dkv: bool):
        self.A.bwd_accumulate(q, k, v, do, prep, dq_acc, dk_acc, dv_acc, causal=causal_flag, scale=scale,
                              first_dq=first_dq, first_dkv=first_dkv)

    def accumulate(self, acc, src, first: bool, out=None):
        self.A.accumulate(acc, src, first=first, out=out)


# ------------------------------------------------------------------ per-rank work
def _check_shards(q, k, v):
    if q.dim() != 5 or k.dim() != 5 or q.shape[0] != 2 or k.shape[0] != 2:
        raise ValueError("shards must be [2, B, H, C, D]")
    if k.shape != v.shape or q.shape[1] != k.shape[1] or q.shape[3:] != k.shape[3:]:
        raise ValueError("q [2,B,Hq,C,D] and k, v [2,B,Hkv,C,D] must agree")


class _Lanes:
    """Two CUDA streams on which the pairs of one ring step that write disjoint
    sums run side by side, so the last, partly filled wave of one pair's
    persistent launch overlaps the start of the other lane's launch.  A step
    runs in rounds; each round forks both lanes from the current stream and
    joins them back into it.  With CPU tensors (the float64 reference ops of
    the tests) the calls simply run in order."""

    def __init__(self, like: torch.Tensor):
        self.streams = [torch.cuda.Stream(like.device), torch.cuda.Stream(like.device)] if like.is_cuda else None

    def run(self, rounds):
        """rounds: [[calls of lane 0, calls of lane 1], ...]"""
        if self.streams is None:
            for rnd in rounds:
                for lane in rnd:
                    for f in lane:
                        f()
            return
        cur = torch.cuda.current_stream(self.streams[0].device)
        for rnd in rounds:
            for st, lane in zip(self.streams, rnd):
                if not lane:
                    continue
                st.wait_stream(cur)
                with torch.cuda.stream(st):
                    for f in lane:
                        f()
            for st, lane in zip(self.streams, rnd):
                if lane:
                    cur.wait_stream(st)


def _last_use(plans) -> dict[int, tuple[int, int]]:
    last = {}
    for s, (_, pairs) in enumerate(plans):
        for i, (qs, _, _) in enumerate(pairs):
            last[qs] = (s, i)
    if set(last) != {0, 1}:
        raise RuntimeError("ring plan leaves a query chunk without keys")
    return last


class _FwdRank:
    """One rank's forward: running (O, LSE) of its two query chunks."""

    def __init__(self, ops, rank, world, q, causal, scale):
        self.ops, self.q, self.scale = ops, q, scale
        self.plans = ring_plans(rank, world, causal)
        self.last = _last_use(self.plans)
        self.o_acc = ops.empty_acc(q.shape, q)
        self.lse = ops.empty_acc(q.shape[:-1], q)
        self.out = torch.empty_like(q)
        self.started = [False, False]
        self.lanes = _Lanes(q)

    def step(self, s, k_cur, v_cur):
        # the pairs of query chunk qs fold into its own running result: lane qs
        lanes = [[], []]
        for i, (qs, ks, cflag) in enumerate(self.plans[s][1]):
            lanes[qs].append(functools.partial(
                self.ops.fwd_merge, self.q[qs], k_cur[ks], v_cur[ks], cflag, self.scale, self.o_acc[qs],
                self.lse[qs], first=not self.started[qs], out=self.out[qs] if self.last[qs] == (s, i) else None))
            self.started[qs] = True
        self.lanes.run([lanes])


class _BwdRank:
    """One rank's backward: row statistics once per query chunk, local fp32
    dQ sums, pair gradients added straight into the travelling dK/dV sums."""

    def __init__(self, ops, rank, world, q, o, do, lse, causal, scale):
        self.ops, self.q, self.do, self.scale = ops, q, do, scale
        # fa_bwd_stats reads LSE one element at a time (4-byte alignment)
        self.prep = [ops.bwd_prepare(o[i], do[i], lse[i], scale) for i in (0, 1)]
        self.plans = ring_plans(rank, world, causal)
        self.last = _last_use(self.plans)
        self.dq_acc = ops.empty_acc(q.shape, q)
        self.dq = torch.empty_like(q)
        self.started = [False, False]
        self.lanes = _Lanes(q)

    def step(self, s, k_cur, v_cur, dk_acc, dv_acc):
        """Step s's pairs: dQ into the local sums, dK/dV into the sums of the
        shard this rank holds (fresh at step 0, when the shard is its own).
        Pair (qs, ks) writes the sums of query chunk qs and key chunk ks, so
        the pairs run in two rounds, (0,0) beside (1,1), then (0,1) beside
        (1,0): lane qs, and no two pairs of a round share a sum.  The first /
        last flags follow that execution order."""
        pairs = self.plans[s][1]
        order = [e for r in (0, 1) for e in enumerate(pairs) if (e[1][0] + e[1][1]) % 2 == r]
        final = {qs: max(pos for pos, (_, (q2, _, _)) in enumerate(order) if q2 == qs)
                 for qs in (0, 1) if self.last[qs][0] == s}
        rounds = [[[], []], [[], []]]
        touched = [False, False]
        for pos, (i, (qs, ks, cflag)) in enumerate(order):
            lane = rounds[(qs + ks) % 2][qs]
            lane.append(functools.partial(
                self.ops.bwd_accumulate, self.q[qs], k_cur[ks], v_cur[ks], self.do[qs], self.prep[qs], cflag,
                self.scale, self.dq_acc[qs], dk_acc[ks], dv_acc[ks], first_dq=not self.started[qs],
                first_dkv=s == 0 and not touched[ks]))
            self.started[qs] = True
            touched[ks] = True
            if final.get(qs) == pos:
                lane.append(functools.partial(self.ops.accumulate, self.dq_acc[qs], None, first=False,
                                              out=self.dq[qs]))
        self.lanes.run(rounds)
        if s == 0:
            for ks in (0, 1):
                if not touched[ks]:
                    self.ops.accumulate(dk_acc[ks], None, first=True)
                    self.ops.accumulate(dv_acc[ks], None, first=True)


def _default_scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


# ------------------------------------------------------------------ all ranks in one process
def virtual_ring_fwd(q_shards, k_shards, v_shards, causal: bool = True, scale: float | None = None, ops=None):
    """The ring forward of len(q_shards) ranks run in one process (one device),
    shard by shard in the ring's own order: the same pairs, merges and
    arithmetic as ring_attention_fwd, with the exchange replaced by indexing.
    Returns [(o shard, lse shard)] per rank."""
    ops = KernelOps() if ops is None else ops
    R = len(q_shards)
    for r in range(R):
        _check_shards(q_shards[r], k_shards[r], v_shards[r])
    scale = _default_scale(q_shards[0], scale)
    ranks = [_FwdRank(ops, r, R, q_shards[r], causal, scale) for r in range(R)]
    for s in range(R):
        for r in range(R):
            src = (r - s) % R
            ranks[r].step(s, k_shards[src], v_shards[src])
    return [(rk.out, rk.lse) for rk in ranks]


def virtual_ring_bwd(q_shards, k_shards, v_shards, o_shards, do_shards, lse_shards, causal: bool = True,
                     scale: float | None = None, ops=None):
    """The ring backward of len(q_shards) ranks in one process; the dK/dV sums
    of shard `src` receive their terms in the same order as on the ring
    (rank src at step 0, rank src+1 at step 1, ...).  Returns [(dq, dk, dv)]."""
    ops = KernelOps() if ops is None else ops
    R = len(q_shards)
    scale = _default_scale(q_shards[0], scale)
    ranks = [_BwdRank(ops, r, R, q_shards[r], o_shards[r], do_shards[r], lse_shards[r], causal, scale)
             for r in range(R)]
    dk_acc = [ops.empty_acc(k.shape, k) for k in k_shards]
    dv_acc = [ops.empty_acc(v.shape, v) for v in v_shards]
    for s in range(R):
        for r in range(R):
            src = (r - s) % R
            ranks[r].step(s, k_shards[src], v_shards[src], dk_acc[src], dv_acc[src])
    out = []
    for r in range(R):
        dk, dv = torch.empty_like(k_shards[r]), torch.empty_like(v_shards[r])
        ops.accumulate(dk_acc[r], None, first=False, out=dk)
        ops.accumulate(dv_acc[r], None, first=False, out=dv)
        out.append((ranks[r].dq, dk, dv))
    return out


# ------------------------------------------------------------------ the ring over torch.distributed
class _RingComm:
    """Send to rank r+1 and receive from rank r-1 of `group` (batched P2P)."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        to_global = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
        self.next = to_global((self.rank + 1) % self.world)
        self.prev = to_global((self.rank - 1) % self.world)

    def shift(self, tensors, into):
        """Post the transfer; returns the works to wait on (send and receive)."""
        p2p = []
        for t, buf in zip(tensors, into):
            p2p.append(dist.P2POp(dist.isend, t, self.next, self.group))
            p2p.append(dist.P2POp(dist.irecv, buf, self.prev, self.group))
        return dist.batch_isend_irecv(p2p)


def _wait(works):
    for w in works:
        w.wait()


def ring_attention_fwd(q, k, v, causal: bool = True, scale: float | None = None, group=None, ops=None):
    """This rank's part of the attention of a zigzag-sharded sequence.

    q [2, B, Hq, C, D], k, v [2, B, Hkv, C, D]: this rank's shards
    (shard_sequence).  Every rank of `group` calls this with its own shards.
    Returns (o [2, B, Hq, C, D], lse [2, B, Hq, C]) of this rank's queries
    over the whole sequence."""
    ops = KernelOps() if ops is None else ops
    _check_shards(q, k, v)
    comm = _RingComm(group)
    R = comm.world
    scale = _default_scale(q, scale)
    me = _FwdRank(ops, comm.rank, R, q, causal, scale)
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2 if R > 2 else min(R - 1, 1))]
    cur = (k, v)
    for s in range(R):
        works = comm.shift(cur, bufs[s % 2]) if s + 1 < R else None
        me.step(s, *cur)
        if works is not None:
            _wait(works)
            cur = bufs[s % 2]
    return me.out, me.lse


def ring_attention_bwd(q, k, v, o, do, lse, causal: bool = True, scale: float | None = None, group=None,
                       ops=None):
    """Gradients of this rank's shards: (dq [2,B,Hq,C,D], dk, dv [2,B,Hkv,C,D]).
    o and lse are this rank's outputs of ring_attention_fwd (the full rows'
    statistics); do is the incoming gradient of o."""
    ops = KernelOps() if ops is None else ops
    _check_shards(q, k, v)
    comm = _RingComm(group)
    R = comm.world
    scale = _default_scale(q, scale)
    me = _BwdRank(ops, comm.rank, R, q, o, do, lse, causal, scale)
    n_kv = 2 if R > 2 else min(R - 1, 1)
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(n_kv)]
    acc = [(ops.empty_acc(k.shape, k), ops.empty_acc(v.shape, v)) for _ in range(2 if R > 1 else 1)]
    cur = (k, v)
    acc_cur = acc[0]
    acc_works = None
    for s in range(R):
        kv_works = comm.shift(cur, kv_bufs[s % 2]) if s + 1 < R else None
        if acc_works is not None:
            _wait(acc_works)
            acc_cur = acc[s % 2]
        me.step(s, *cur, *acc_cur)
        if R > 1:
            # the sums move on every step, the last hop bringing them home
            acc_works = comm.shift(acc_cur, acc[(s + 1) % 2])
        if kv_works is not None:
            _wait(kv_works)
            cur = kv_bufs[s % 2]
    if acc_works is not None:
        _wait(acc_works)
        acc_cur = acc[R % 2]
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    ops.accumulate(acc_cur[0], None, first=False, out=dk)
    ops.accumulate(acc_cur[1], None, first=False, out=dv)
    return me.dq, dk, dv
