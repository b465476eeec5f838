"""The fused steps of sequence-sharded attention against the fp64 oracle.

fa_fwd_merge folds one key block's attention into a running fp32 result in
the forward kernel's epilogue; fa_bwd_stats + fa_bwd_accumulate form a query
block's row statistics once and add each key block's gradient terms into fp32
sums in the backward kernels' epilogues.  Here a query block of N rows meets
two key blocks of N keys each (the first "below the diagonal": unmasked, the
second "on it": causal), exactly the pairs a context-parallel rank computes,
and the merged / summed results are compared with the oracle's block
functions joined by its log-sum-exp merge (oracle.attention_forward_block,
merge_partials, attention_backward_block), at the parity tolerances.  The
backward steps run in both backward modes: the fused kernel (default for
D = 128; dQ reduced straight into the fp32 sum) and the separate passes.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, G_TOL = 2e-2, 1e-3, 2e-2


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * math.sqrt(b.size)))


def _f64(t):
    return t.float().cpu().double().numpy()


@pytest.mark.parametrize("mode", ["auto", "deterministic"])
@pytest.mark.parametrize("B,Hq,Hkv,N,D", [(1, 4, 2, 300, 128), (2, 2, 2, 256, 64), (1, 8, 1, 1000, 128)])
def test_fused_pair_steps_match_oracle(B, Hq, Hkv, N, D, mode):
    dev = _gpu()
    with A.bwd_mode(mode):
        _pair_steps(dev, B, Hq, Hkv, N, D)


def _pair_steps(dev, B, Hq, Hkv, N, D):
    g = torch.Generator().manual_seed(4000 + N + D)
    q, do = (torch.randn(B, Hq, N, D, generator=g).to(torch.bfloat16) for _ in range(2))
    k0, v0, k1, v1 = (torch.randn(B, Hkv, N, D, generator=g).to(torch.bfloat16) for _ in range(4))
    sc = 1.0 / math.sqrt(D)
    # oracle: the query block sits at offset N, key block 0 at 0 (unmasked), key block 1 at N (diagonal)
    o0, l0 = oracle.attention_forward_block(q, k0, v0, sc, True, N, 0)
    o1, l1 = oracle.attention_forward_block(q, k1, v1, sc, True, N, N)
    o_ref, lse_ref = oracle.merge_partials([o0, o1], [l0, l1])

    qd, dod, k0d, v0d, k1d, v1d = (x.to(dev) for x in (q, do, k0, v0, k1, v1))
    o_acc = torch.empty(B, Hq, N, D, device=dev, dtype=torch.float32)
    lse_acc = torch.empty(B, Hq, N, device=dev, dtype=torch.float32)
    out = torch.empty(B, Hq, N, D, device=dev, dtype=torch.bfloat16)
    A.fwd_merge(qd, k0d, v0d, o_acc, lse_acc, causal=False, scale=sc, first=True)
    A.fwd_merge(qd, k1d, v1d, o_acc, lse_acc, causal=True, scale=sc, first=False, out=out)
    assert A.device_status(dev) == A.FA_OK
    assert np.abs(_f64(o_acc) - o_ref).max() <= O_TOL
    assert np.abs(_f64(out) - o_ref).max() <= O_TOL
    assert np.abs(_f64(lse_acc) - lse_ref).max() <= LSE_TOL

    # backward of the same pairs: statistics of the query block once, two accumulating calls
    dq0, dk0, dv0 = oracle.attention_backward_block(q, k0, v0, o_ref, do, lse_ref, sc, True, N, 0)
    dq1, dk1, dv1 = oracle.attention_backward_block(q, k1, v1, o_ref, do, lse_ref, sc, True, N, N)
    ws = A.bwd_stats(out, dod, lse_acc, scale=sc)
    dq_acc = torch.full((B, Hq, N, D), float("nan"), device=dev)      # overwritten by the first call
    dk_acc = [torch.full((B, Hkv, N, D), float("nan"), device=dev) for _ in range(2)]
    dv_acc = [torch.full((B, Hkv, N, D), float("nan"), device=dev) for _ in range(2)]
    A.bwd_accumulate(qd, k0d, v0d, dod, ws, dq_acc, dk_acc[0], dv_acc[0], causal=False, scale=sc,
                     first_dq=True, first_dkv=True)
    A.bwd_accumulate(qd, k1d, v1d, dod, ws, dq_acc, dk_acc[1], dv_acc[1], causal=True, scale=sc,
                     first_dq=False, first_dkv=True)
    # adding (not first) into existing sums: a second pass over block 0 doubles its terms
    A.bwd_accumulate(qd, k0d, v0d, dod, ws, dq_acc, dk_acc[0], dv_acc[0], causal=False, scale=sc,
                     first_dq=False, first_dkv=False)
    assert A.device_status(dev) == A.FA_OK
    for name, got, ref in (("dq", dq_acc, 2 * dq0 + dq1), ("dk0", dk_acc[0], 2 * dk0), ("dv0", dv_acc[0], 2 * dv0),
                           ("dk1", dk_acc[1], dk1), ("dv1", dv_acc[1], dv1)):
        e = rel_fro(_f64(got), ref)
        assert e <= G_TOL, f"{name} rel err {e}"
