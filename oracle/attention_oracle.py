"""fp64 CPU oracle for exact (tiled) scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library and imports nothing from it; the product path never
calls it.

Everything here is computed in float64 from the exact bf16 input values.  The
functions are the plain definitions, written so that they can be checked
against the pages by eye:

* Standard attention (FlashAttention V2 deep dive, section "Attention反向传播的
  「内存泄漏」难题", the standard-forward listing; Ascend ops-transformer
  article, section 一 "标准注意力"):  S = Q K^T * scale, P = softmax(S) row-wise,
  O = P V.  The per-row log-sum-exp  lse_i = log sum_j exp(s_ij)  is the
  statistic the forward hands to the backward (deep dive, section 改进3,
  "log-sum-exp 的计算顺序").
* Backward by recomputation (deep dive, section 改进1 "IO感知的算子调度"):
  P is recomputed from the saved statistic instead of being stored.  The
  gradient of the softmax is the closed form  dS = P o (dP - D),
  D_i = sum_j P_ij dP_ij.  The listing on that page multiplies dP by
  (P - P^2), which is only the diagonal of the softmax Jacobian; the closed
  form is used instead (the listing's rule is kept as a negative test).
* The blocked variant (FlashAttention glossary, sections 2.1 "分块计算", 2.2
  "在线Softmax", 2.3 "完整算法流程"; Ascend article, section 三 "增量 Softmax"):
  Q is cut into row blocks, K/V into column blocks, and a running max m and
  running sum l per row are updated block by block with the final O / l
  correction.  The glossary's listing leaves the inner loop over j implicit,
  takes the block max over all rows at once, and rescales O by a factor that
  is always 1; this variant follows the per-row update the prose describes.

Conventions: q, do are [B, Hq, N, D]; k, v are [B, Hkv, N, D]; query head h
reads K/V head h // (Hq // Hkv) (contiguous groups).  Causal means key j is
visible to query i iff j <= i (for Nq new queries over an Nk-long K/V
history, attention_forward_kv: iff j <= Nk - Nq + i).  lse is the natural log
of the scaled logits.
Parity status: every function here is pinned, by tests/test_oracle_pins.py
(closed forms, invariants, hand-worked golden values, brute force, central
finite differences and a torch autograd cross-check) and, for the
sequence-sharded pieces at the end, tests/test_oracle_sequence_shards.py
(a hand-worked merge, scalar brute force, key and query partitions against
the full-sequence functions above, and a planted mistake).
"""
from __future__ import annotations

import numpy as np

_ROW_CHUNK = 256


def kv_head_of(hq: int, Hq: int, Hkv: int) -> int:
    """GQA head map: contiguous groups of Hq/Hkv query heads share a K/V head."""
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return hq // (Hq // Hkv)


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (possibly bf16)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def scores(q_rows: np.ndarray, k: np.ndarray, scale: float, rows: np.ndarray, causal: bool) -> np.ndarray:
    """s_ij = scale * q_i . k_j for the given query rows; -inf where j > i (causal)."""
    s = scale * (q_rows @ k.T)
    if causal:
        cols = np.arange(k.shape[0])
        s = np.where(cols[None, :] > rows[:, None], -np.inf, s)
    return s


def row_lse(s: np.ndarray) -> np.ndarray:
    """lse_i = log sum_j exp(s_ij), evaluated as m_i + log sum_j exp(s_ij - m_i)."""
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


def probs(s: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """p_ij = exp(s_ij - lse_i)  (row-wise softmax of the scaled logits)."""
    return np.exp(s - lse[:, None])


def _head_forward(qh, kh, vh, scale, causal, rows=None):
    N = kh.shape[0]
    rows = np.arange(qh.shape[0]) if rows is None else np.asarray(rows)
    o = np.empty((len(rows), vh.shape[1]))
    lse = np.empty(len(rows))
    for c0 in range(0, len(rows), _ROW_CHUNK):
        r = rows[c0:c0 + _ROW_CHUNK]
        s = scores(qh[r], kh, scale, r, causal)
        l = row_lse(s)
        p = probs(s, l)
        o[c0:c0 + len(r)] = p @ vh
        lse[c0:c0 + len(r)] = l
    assert N == kh.shape[0]
    return o, lse


def attention_forward(q, k, v, scale: float, causal: bool):
    """Naive attention, every (b, h): returns (O [B,Hq,N,D], LSE [B,Hq,N]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            o[b, h], lse[b, h] = _head_forward(q[b, h], k[b, g], v[b, g], scale, causal)
    return o, lse


def attention_forward_kv(q, k, v, scale: float, causal: bool):
    """Attention of Nq new queries over an Nk-long K/V history (Nq <= Nk).

    This is the incremental computation with a reused KV cache that the
    Ascend ops-transformer article lists among FlashAttention's suitable cases
    (section 七, multi-turn dialogue).  The pages fix no mask convention for
    it; the plainest reading is used: the new queries are the last Nq
    positions of the sequence, so query i stands at position Nk - Nq + i and,
    with causal masking, sees keys j <= Nk - Nq + i.  With Nq == Nk this is
    attention_forward.  q [B, Hq, Nq, D]; k, v [B, Hkv, Nk, D].  Returns
    (O [B, Hq, Nq, D], LSE [B, Hq, Nq]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    if Nq > Nk:
        raise ValueError("need Nq <= Nk")
    pos = np.arange(Nq) + (Nk - Nq)  # absolute positions of the queries
    o = np.empty_like(q)
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for c0 in range(0, Nq, _ROW_CHUNK):
                sl = slice(c0, min(Nq, c0 + _ROW_CHUNK))
                s = scores(q[b, h, sl], k[b, g], scale, pos[sl], causal)
                l = row_lse(s)
                o[b, h, sl] = probs(s, l) @ v[b, g]
                lse[b, h, sl] = l
    return o, lse


def attention_forward_rows(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """O and LSE of the listed query rows of head (b, h) only (same definition)."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = kv_head_of(h, Hq, Hkv)
    return _head_forward(_f64(q[b, h]), _f64(k[b, g]), _f64(v[b, g]), scale, causal, rows)


def _head_backward(qh, kh, vh, doh, scale, causal, dk_acc, dv_acc, rows=None):
    """Closed-form gradients of L = <O, dO> for one query head.

    dV_j += sum_i p_ij dO_i;  dP_ij = dO_i . v_j;  D_i = sum_j p_ij dP_ij;
    dS_ij = p_ij (dP_ij - D_i);  dQ_i = scale sum_j dS_ij k_j;
    dK_j += scale sum_i dS_ij q_i.
    With `rows` given, only those query rows contribute (their dQ rows are
    returned, in order, and their terms are added to dK/dV); by default all.
    """
    rows = np.arange(qh.shape[0]) if rows is None else np.asarray(rows)
    dq = np.empty((len(rows), qh.shape[1]))
    for c0 in range(0, len(rows), _ROW_CHUNK):
        r = rows[c0:c0 + _ROW_CHUNK]
        s = scores(qh[r], kh, scale, r, causal)
        p = probs(s, row_lse(s))
        dp = doh[r] @ vh.T
        Di = (p * dp).sum(axis=1)
        ds = p * (dp - Di[:, None])
        dq[c0:c0 + len(r)] = scale * (ds @ kh)
        dk_acc += scale * (ds.T @ qh[r])
        dv_acc += p.T @ doh[r]
    return dq


def attention_backward(q, k, v, do, scale: float, causal: bool):
    """Gradients (dQ, dK, dV) of L = <Attention(Q,K,V), dO>, fp64.

    GQA: dK/dV of a K/V head are summed over the query heads of its group.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            dq[b, h] = _head_backward(q[b, h], k[b, g], v[b, g], do[b, h], scale, causal, dk[b, g], dv[b, g])
    return dq, dk, dv


def attention_rows_fwd_bwd(q, k, v, do, scale: float, causal: bool, b: int, h: int, rows):
    """Forward and backward terms of the listed query rows of head (b, h):
    (o_rows, lse_rows, dq_rows, dk_part, dv_part), where dk_part/dv_part are
    the contributions of those rows to dK/dV of the head's K/V head.  Summing
    the parts over a partition of the rows gives the full dK/dV."""
    Hq, Hkv = q.shape[1], k.shape[1]
    g = kv_head_of(h, Hq, Hkv)
    qh, kh, vh, doh = _f64(q[b, h]), _f64(k[b, g]), _f64(v[b, g]), _f64(do[b, h])
    o_r, lse_r = _head_forward(qh, kh, vh, scale, causal, rows)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    dq_r = _head_backward(qh, kh, vh, doh, scale, causal, dk, dv, rows)
    return o_r, lse_r, dq_r, dk, dv


def head_row_stats(qh, kh, vh, doh, scale: float, causal: bool):
    """Per-row (lse_i, D_i) of one query head, every row, with D_i = sum_j p_ij dP_ij."""
    N = qh.shape[0]
    lse = np.empty(N)
    Dv = np.empty(N)
    for c0 in range(0, N, _ROW_CHUNK):
        r = np.arange(c0, min(N, c0 + _ROW_CHUNK))
        kcols = (r[-1] + 1) if causal else kh.shape[0]  # columns past the last row are masked anyway
        s = scores(qh[r], kh[:kcols], scale, r, causal)
        l = row_lse(s)
        p = probs(s, l)
        dp = doh[r] @ vh[:kcols].T
        lse[r] = l
        Dv[r] = (p * dp).sum(axis=1)
    return lse, Dv


def attention_backward_sampled(q, k, v, do, scale: float, causal: bool, b: int, hkv: int, q_rows, kv_rows):
    """Sampled gradients for K/V head (b, hkv) and its query-head group.

    Returns (dq [G, len(q_rows), D], dk [len(kv_rows), D], dv [len(kv_rows), D]),
    where G = Hq/Hkv query heads of the group in order.  Column j of the
    gradient needs p_ij and D_i for every row i, so the full per-row
    statistics of each head are computed first (head_row_stats).
    """
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    kh, vh = _f64(k[b, hkv]), _f64(v[b, hkv])
    q_rows = np.asarray(q_rows)
    kv_rows = np.asarray(kv_rows)
    N = kh.shape[0]
    dq = np.empty((G, len(q_rows), kh.shape[1]))
    dk = np.zeros((len(kv_rows), kh.shape[1]))
    dv = np.zeros((len(kv_rows), kh.shape[1]))
    for gi in range(G):
        h = hkv * G + gi
        qh, doh = _f64(q[b, h]), _f64(do[b, h])
        lse, Dv = head_row_stats(qh, kh, vh, doh, scale, causal)
        # dQ rows: dQ_i = scale * sum_j p_ij (dP_ij - D_i) k_j
        s = scores(qh[q_rows], kh, scale, q_rows, causal)
        p = probs(s, lse[q_rows])
        dp = doh[q_rows] @ vh.T
        dq[gi] = scale * ((p * (dp - Dv[q_rows][:, None])) @ kh)
        # dK/dV columns: need every row i (all rows i >= j when causal)
        allr = np.arange(N)
        sc = scale * (qh @ kh[kv_rows].T)  # [N, J]
        if causal:
            sc = np.where(kv_rows[None, :] > allr[:, None], -np.inf, sc)
        pc = np.exp(sc - lse[:, None])
        dpc = doh @ vh[kv_rows].T
        dsc = pc * (dpc - Dv[:, None])
        dk += scale * (dsc.T @ qh)
        dv += pc.T @ doh
    return dq, dk, dv


def attention_forward_blocked(q, k, v, scale: float, causal: bool, block_r: int = 64, block_c: int = 64):
    """Tiled forward with the online (incremental) softmax, fp64.

    For each row block Q_i and each column block K_j, V_j:
      S_ij = scale Q_i K_j^T (masked);  m_new = max(m, rowmax S_ij);
      P~ = exp(S_ij - m_new);  l = exp(m - m_new) l + rowsum P~;
      O = exp(m - m_new) O + P~ V_j;  m = m_new.
    Finally O = O / l and lse = m + log l.  Block sizes need not divide N.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            kh, vh = k[b, g], v[b, g]
            for i0 in range(0, N, block_r):
                rows = np.arange(i0, min(N, i0 + block_r))
                qi = q[b, h, rows]
                m = np.full(len(rows), -np.inf)
                l = np.zeros(len(rows))
                acc = np.zeros((len(rows), D))
                for j0 in range(0, N, block_c):
                    cols = np.arange(j0, min(N, j0 + block_c))
                    if causal and cols[0] > rows[-1]:
                        break  # block entirely above the diagonal
                    s = scale * (qi @ kh[cols].T)
                    if causal:
                        s = np.where(cols[None, :] > rows[:, None], -np.inf, s)
                    m_new = np.maximum(m, s.max(axis=1))
                    pt = np.exp(s - m_new[:, None])
                    alpha = np.exp(m - m_new)
                    l = alpha * l + pt.sum(axis=1)
                    acc = alpha[:, None] * acc + pt @ vh[cols]
                    m = m_new
                o[b, h, rows] = acc / l[:, None]
                lse[b, h, rows] = m + np.log(l)
    return o, lse


# ---------------------------------------------------------------------------
# Sequence-sharded attention (FlashAttention glossary, section 3.2 "FlashAttention
# v2改进", item 2 "序列并行"): the sequence is split across devices and each
# device works on its part.  The page says the per-device attention results
# are summed (AllReduce); a plain sum of the per-shard outputs is not the
# attention of the whole sequence.  What is exact is the log-sum-exp merge
# below: a shard's result over a block of keys is the softmax restricted to
# those keys, and re-weighting each by the share of the row's total exp-mass
# that falls in its block gives the full softmax.  The functions here are that
# definition written out for one key block at a time; positions are absolute
# (q_off, k_off), so causal masking compares the rows' and keys' places in the
# whole sequence.


def _block_mask(n_q: int, n_k: int, q_off: int, k_off: int, causal: bool) -> np.ndarray:
    """visible[i, j]: key k_off + j may be seen by query q_off + i."""
    if not causal:
        return np.ones((n_q, n_k), dtype=bool)
    return (np.arange(n_k)[None, :] + k_off) <= (np.arange(n_q)[:, None] + q_off)


def attention_forward_block(q, k, v, scale: float, causal: bool, q_off: int = 0, k_off: int = 0):
    """Attention of the queries q (absolute positions q_off ...) over ONE block
    of keys k, v (positions k_off ...), normalised over that block only.

    Returns (O_part [B,Hq,Nq,D], LSE_part [B,Hq,Nq]) in fp64 with
    LSE_part_i = log sum_{j in block, visible} exp(s_ij) and
    O_part_i = sum_j exp(s_ij - LSE_part_i) v_j.  A row that sees no key of
    the block gets O_part = 0 and LSE_part = -inf (it carries no mass)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    vis = _block_mask(Nq, Nk, q_off, k_off, causal)
    o = np.zeros_like(q)
    lse = np.full((B, Hq, Nq), -np.inf)
    seen = vis.any(axis=1)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            for c0 in range(0, Nq, _ROW_CHUNK):
                sl = slice(c0, min(Nq, c0 + _ROW_CHUNK))
                rows = np.nonzero(seen[sl])[0] + c0
                if len(rows) == 0:
                    continue
                s = scale * (q[b, h, rows] @ k[b, g].T)
                s = np.where(vis[rows], s, -np.inf)
                l = row_lse(s)
                o[b, h, rows] = probs(s, l) @ v[b, g]
                lse[b, h, rows] = l
    return o, lse


def merge_partials(o_parts, lse_parts):
    """Combine the partial results of disjoint key blocks into the result over
    their union:  LSE = log sum_r exp(LSE_r),  O = sum_r exp(LSE_r - LSE) O_r.

    o_parts: sequence of [..., D] arrays; lse_parts: matching [...] arrays.
    Rows whose every part is -inf stay O = 0, LSE = -inf."""
    lse_stack = np.stack([_f64(x) for x in lse_parts])
    o_stack = np.stack([_f64(x) for x in o_parts])
    m = lse_stack.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w_raw = np.exp(lse_stack - m_safe[None])          # 0 for -inf parts
    total = w_raw.sum(axis=0)
    lse = np.where(total > 0, m_safe + np.log(np.where(total > 0, total, 1.0)), -np.inf)
    w = np.where(total[None] > 0, w_raw / np.where(total > 0, total, 1.0)[None], 0.0)
    o = (w[..., None] * o_stack).sum(axis=0)
    return o, lse


def attention_backward_block(q, k, v, o, do, lse, scale: float, causal: bool, q_off: int = 0, k_off: int = 0):
    """Gradient terms of L = <O, dO> that involve ONE block of keys, given the
    whole rows' statistics: o (the full attention output) and lse (the full
    log-sum-exp), as the recomputation of the deep dive's section 改进1 uses
    them.  With p_ij = exp(s_ij - lse_i) over the block's visible keys:
        dV_j = sum_i p_ij dO_i,   dP_ij = dO_i . v_j,   D_i = dO_i . o_i,
        dS_ij = p_ij (dP_ij - D_i),
        dQ_i^(block) = scale sum_{j in block} dS_ij k_j,   dK_j = scale sum_i dS_ij q_i.
    D_i = dO_i . o_i equals sum over ALL keys of p_ij dP_ij because
    o_i = sum_j p_ij v_j.  Summing dQ^(block) over a partition of the keys gives
    dQ; dK, dV of a key come from its own block alone (summed over the query
    blocks and over a GQA group's query heads).
    Returns (dQ_part [B,Hq,Nq,D], dK [B,Hkv,Nk,D], dV [B,Hkv,Nk,D]) in fp64."""
    q, k, v, o, do, lse = _f64(q), _f64(k), _f64(v), _f64(o), _f64(do), _f64(lse)
    B, Hq, Nq, D = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    vis = _block_mask(Nq, Nk, q_off, k_off, causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            kh, vh = k[b, g], v[b, g]
            for c0 in range(0, Nq, _ROW_CHUNK):
                r = np.arange(c0, min(Nq, c0 + _ROW_CHUNK))
                s = np.where(vis[r], scale * (q[b, h, r] @ kh.T), -np.inf)
                p = np.exp(s - lse[b, h, r][:, None])
                dp = do[b, h, r] @ vh.T
                Di = (do[b, h, r] * o[b, h, r]).sum(axis=1)
                ds = p * (dp - Di[:, None])
                dq[b, h, r] = scale * (ds @ kh)
                dk[b, g] += scale * (ds.T @ q[b, h, r])
                dv[b, g] += p.T @ do[b, h, r]
    return dq, dk, dv
