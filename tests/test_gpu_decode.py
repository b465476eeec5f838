"""GPU parity of fa_decode (Nq new queries over an Nk-long K/V history,
split over the key axis) against the fp64 oracle's attention_forward_kv.

Inputs are bf16 and the kernel rounds P to bf16 for the P V product, as the
square forward does, so the forward tolerances apply:
  O max abs <= 2e-2, LSE max abs <= 1e-3.
Shapes cover one and several key ranges, partial last key tiles, GQA groups
whose rows span several 16-row blocks, Nq == Nk, both masks and D = 64, 128.
"""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import KV_WORKLOADS, KvWorkload, make_kv_inputs

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-3


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


SMALL = [
    # B, Hq, Hkv, Nq, Nk, D, causal
    (1, 2, 2, 1, 1, 128, True),
    (1, 2, 2, 1, 200, 128, True),
    (2, 8, 2, 1, 1000, 128, True),
    (1, 8, 1, 3, 777, 64, True),      # 24 rows per K/V head: two row blocks
    (1, 4, 4, 16, 100, 128, True),
    (1, 2, 2, 5, 5, 128, True),       # Nq == Nk: the square causal case
    (1, 16, 2, 2, 4096, 128, False),
    (1, 2, 1, 17, 300, 64, True),
    (3, 4, 2, 4, 9000, 128, True),    # many key ranges
    (1, 64, 8, 1, 129, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,D,causal", SMALL)
def test_decode_small(B, Hq, Hkv, Nq, Nk, D, causal):
    dev = _gpu()
    wl = KvWorkload("dec", B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, D=D, causal=causal, seed=3000 + Nk + Nq)
    q, k, v = make_kv_inputs(wl)
    o, lse = A.decode(q.to(dev), k.to(dev), v.to(dev), causal=causal)
    assert A.device_status(dev) == A.FA_OK, f"sites {A.timeout_sites():#x}"
    o_ref, lse_ref = oracle.attention_forward_kv(q, k, v, wl.softmax_scale, causal)
    eo = np.abs(o.float().cpu().double().numpy() - o_ref).max()
    el = np.abs(lse.double().cpu().numpy() - lse_ref).max()
    assert eo <= O_TOL, f"O max abs err {eo}"
    assert el <= LSE_TOL, f"LSE max abs err {el}"


def test_decode_matches_last_rows_of_square_kernel():
    """The suffix identity on the GPU: decoding the last Nq queries equals the
    last Nq rows of the square causal forward kernel (two independent
    kernels; bf16 outputs compared at the parity tolerance)."""
    dev = _gpu()
    wl = KvWorkload("suffix", B=1, Hq=8, Hkv=2, Nq=1000, Nk=1000, D=128, causal=True, seed=41)
    q, k, v = (x.to(dev) for x in make_kv_inputs(wl))
    o_sq, lse_sq = A.fwd(q, k, v, causal=True)
    for nq in (1, 7, 64):
        o, lse = A.decode(q[:, :, -nq:].contiguous(), k, v, causal=True)
        assert (o.float() - o_sq[:, :, -nq:].float()).abs().max().item() <= O_TOL
        assert (lse - lse_sq[:, :, -nq:]).abs().max().item() <= LSE_TOL


@pytest.mark.timeout(900)
def test_decode_workload_full_size():
    """The bench configuration (B=8, 64 query over 8 K/V heads, Nk=32768),
    launched in full; every query row of three (batch, K/V head) groups
    checked against the oracle, the rest for finiteness."""
    dev = _gpu()
    wl = KV_WORKLOADS["decode70b"]
    q, k, v = make_kv_inputs(wl)
    o, lse = A.decode(q.to(dev), k.to(dev), v.to(dev), causal=wl.causal)
    assert A.device_status(dev) == A.FA_OK
    o = o.float().cpu().double().numpy()
    lse = lse.double().cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    G = wl.Hq // wl.Hkv
    for b, hk in ((0, 0), (3, 5), (7, 7)):
        hs = slice(hk * G, (hk + 1) * G)
        o_ref, lse_ref = oracle.attention_forward_kv(q[b:b + 1, hs], k[b:b + 1, hk:hk + 1], v[b:b + 1, hk:hk + 1],
                                                     wl.softmax_scale, wl.causal)
        assert np.abs(o[b, hs] - o_ref[0]).max() <= O_TOL
        assert np.abs(lse[b, hs] - lse_ref[0]).max() <= LSE_TOL


def test_decode_repeat_calls_identical():
    """No reductions with varying order: repeated calls are bitwise equal."""
    dev = _gpu()
    wl = KvWorkload("rep", B=2, Hq=8, Hkv=2, Nq=2, Nk=5000, D=128, causal=True, seed=9)
    q, k, v = (x.to(dev) for x in make_kv_inputs(wl))
    a = A.decode(q, k, v)
    b = A.decode(q, k, v)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
