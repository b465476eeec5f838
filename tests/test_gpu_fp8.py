"""GPU parity of the FP8 (e4m3) forward against the fp64 oracle.

The oracle is the plain attention definition applied to the values the e4m3
tensors stand for (element x descale, widened exactly to fp64); nothing about
FP8 enters its arithmetic.  The kernel differs from that exact result in one
deliberate step: the probabilities P (fp32, <= 2^8 with the kernel's stale
row max) are rounded to e4m3 for the P V product.  Rounding to a 3-bit
mantissa has relative error at most 2^-4 and RMS at most 2^-4 / sqrt(3)
(about 0.036) over a binade; those errors are independent across keys, so the
relative Frobenius error of O is about that RMS whatever the attention
spread.  Tolerances:

  LSE  max abs                      <= 1e-3   (row sums use unrounded fp32 P)
  O    ||O - O_ref||_F / ||O_ref||_F <= 5e-2   (the RMS above, with margin)
  O    max abs                      <= 2^-4 * max|V| + 2^-7
"""

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import WORKLOADS, Workload, make_fp8_inputs

pytestmark = pytest.mark.gpu

LSE_TOL, O_REL_TOL = 1e-3, 5e-2


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _dequant(x8, s):
    return x8.to(torch.float64) * s


def _check(o, lse, o_ref, lse_ref, vmax, what):
    el = float(np.abs(lse - lse_ref).max())
    eo = float(np.abs(o - o_ref).max())
    rel = float(np.linalg.norm(o - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert el <= LSE_TOL, f"{what}: LSE max abs err {el}"
    assert rel <= O_REL_TOL, f"{what}: O rel Frobenius err {rel}"
    assert eo <= 2.0 ** -4 * vmax + 2.0 ** -7, f"{what}: O max abs err {eo} (max|V| {vmax})"
    return rel


SMALL = [
    # B, Hq, Hkv, N, causal, sigma_qk
    (1, 2, 2, 128, False, 1.0),
    (1, 2, 2, 128, True, 1.0),
    (2, 3, 3, 17, True, 1.0),
    (1, 4, 2, 300, True, 1.0),
    (1, 2, 2, 1, True, 1.0),
    (1, 2, 2, 1000, False, 1.0),
    (1, 2, 2, 640, True, 3.0),
    (1, 8, 1, 513, True, 1.0),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,sqk", SMALL)
def test_fp8_forward_small(B, Hq, Hkv, N, causal, sqk):
    dev = _gpu()
    wl = Workload("fp8", B=B, Hq=Hq, Hkv=Hkv, N=N, D=128, causal=causal, seed=2000 + N, sigma_qk=sqk)
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(wl)
    sc = wl.softmax_scale
    o, lse = A.fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qs, ks, vs, causal=causal, scale=sc)
    assert A.device_status(dev) == A.FA_OK
    v_deq = _dequant(v8, vs)
    o_ref, lse_ref = oracle.attention_forward(_dequant(q8, qs), _dequant(k8, ks), v_deq, sc, causal)
    _check(o.float().cpu().double().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref,
           float(v_deq.abs().max()), f"{wl}")


@pytest.mark.timeout(900)
@pytest.mark.parametrize("name,heads", [("long", [(0, 0), (1, 31)]), ("llama7b", [(0, 0), (7, 31)]),
                                        ("gqa70b", [(0, 0)])])
def test_fp8_forward_workloads(name, heads):
    """Full-size launch (the configuration bench.py times); all rows of the
    listed (batch, K/V head) groups checked."""
    dev = _gpu()
    wl = WORKLOADS[name]
    q8, k8, v8, qs, ks, vs = make_fp8_inputs(wl)
    sc = wl.softmax_scale
    o, lse = A.fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), qs, ks, vs, causal=wl.causal, scale=sc)
    assert A.device_status(dev) == A.FA_OK
    o = o.float().cpu().double().numpy()
    lse = lse.double().cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    G = wl.Hq // wl.Hkv
    for b, hk in heads:
        hs = slice(hk * G, (hk + 1) * G)
        v_deq = _dequant(v8[b:b + 1, hk:hk + 1], vs)
        o_ref, lse_ref = oracle.attention_forward(_dequant(q8[b:b + 1, hs], qs), _dequant(k8[b:b + 1, hk:hk + 1], ks),
                                                  v_deq, sc, wl.causal)
        _check(o[b, hs], lse[b, hs], o_ref[0], lse_ref[0], float(v_deq.abs().max()), f"{name} b={b} hkv={hk}")


def test_fp8_matches_bf16_kernel_on_exact_values():
    """With power-of-two descales every value the e4m3 tensors stand for is
    also exact in bf16, so both kernels see identical inputs: LSE agrees to
    fp32 accumulation order and O differs only by the e4m3 rounding of P."""
    dev = _gpu()
    wl = Workload("fp8x", B=1, Hq=4, Hkv=4, N=384, D=128, causal=True, seed=77)
    q8, k8, v8, _, _, _ = make_fp8_inputs(wl)
    s2 = 2.0 ** -6
    q, k, v = (_dequant(x, s2).to(torch.bfloat16) for x in (q8, k8, v8))
    assert all(torch.equal(_dequant(x8, s2), x.double()) for x8, x in ((q8, q), (k8, k), (v8, v)))
    o16, lse16 = A.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    o8, lse8 = A.fwd_fp8(q8.to(dev), k8.to(dev), v8.to(dev), s2, s2, s2, causal=True)
    assert A.device_status(dev) == A.FA_OK
    d_lse = (lse16 - lse8).abs().max().item()
    rel = ((o16.float() - o8.float()).norm() / o16.float().norm()).item()
    assert d_lse <= 1e-3, d_lse
    assert rel <= O_REL_TOL, rel
