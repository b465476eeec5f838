"""GPU parity of sequence-sharded (context-parallel) attention.

* fa_lse_merge against the oracle's log-sum-exp merge (fp32 arithmetic:
  1e-5 absolute on O and LSE; the bf16 copy within bf16 rounding), including
  rows with no mass on one or both sides and the `first` form;
* fa_accumulate bit for bit against IEEE fp32 addition done by numpy and the
  round-to-nearest-even bf16 conversion of torch on CPU;
* the ring of R ranks run on one GPU (virtual ranks: the same pairs, kernels,
  merges and accumulations as on R GPUs, the exchange replaced by indexing)
  against the full-sequence oracle at the tolerances of the single-kernel
  path: O max abs <= 2e-2, LSE <= 1e-3, gradients rel Frobenius <= 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200 import context_parallel as cp
from tiled_attention_16_b200.workloads import sample_indices

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, G_TOL = 2e-2, 1e-3, 2e-2


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * math.sqrt(b.size)))


def _f64(t):
    return t.detach().float().cpu().double().numpy()


@pytest.mark.parametrize("D", [64, 128])
def test_lse_merge_kernel(D):
    dev = _gpu()
    g = torch.Generator().manual_seed(40 + D)
    shape = (2, 3, 333)
    o_part = (torch.randn(*shape, D, generator=g) * 2).to(torch.bfloat16)
    o_acc = torch.randn(*shape, D, generator=g, dtype=torch.float32)
    lse_part = torch.randn(*shape, generator=g) * 5
    lse_acc = torch.randn(*shape, generator=g) * 5
    lse_part.view(-1)[::7] = -math.inf      # the part saw no key
    lse_acc.view(-1)[::11] = -math.inf      # nothing merged so far has mass
    lse_part.view(-1)[::77] = -math.inf     # (some rows: neither)
    lse_acc.view(-1)[::77] = -math.inf
    o_ref, lse_ref = oracle.merge_partials([o_acc.double().numpy(), o_part.double().numpy()],
                                           [lse_acc.double().numpy(), lse_part.double().numpy()])
    oa, la = o_acc.to(dev), lse_acc.to(dev)
    out = torch.empty_like(o_part, device=dev)
    A.lse_merge(oa, la, o_part.to(dev), lse_part.to(dev), first=False, out=out)
    assert A.device_status() == A.FA_OK
    la_c = la.cpu().double().numpy()
    assert np.array_equal(np.isneginf(la_c), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    assert np.abs(la_c[fin] - lse_ref[fin]).max() <= 1e-5
    assert np.abs(_f64(oa) - o_ref).max() <= 1e-5
    assert np.abs(_f64(out) - o_ref).max() <= 2.0 ** -8 * np.abs(o_ref).max() + 1e-5
    # first: the running result is set from the part (no-mass rows become 0)
    oa2, la2 = torch.full_like(oa, float("nan")), torch.full_like(la, float("nan"))
    A.lse_merge(oa2, la2, o_part.to(dev), lse_part.to(dev), first=True)
    keep = torch.isfinite(lse_part)[..., None]
    assert torch.equal(oa2.cpu(), torch.where(keep, o_part.float(), torch.zeros(())))
    assert torch.equal(la2.cpu(), lse_part)
    # nothing to merge: no launch, no error
    A.lse_merge(oa[:0], la[:0], o_part.to(dev)[:0], lse_part.to(dev)[:0])


def test_accumulate_kernel_bit_exact():
    dev = _gpu()
    g = torch.Generator().manual_seed(50)
    n = 8 * 12345
    acc = torch.randn(n, generator=g, dtype=torch.float32)
    src = torch.randn(n, generator=g).to(torch.bfloat16)
    want = (acc.numpy() + src.float().numpy()).astype(np.float32)     # IEEE fp32 round-to-nearest adds
    a = acc.to(dev)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    A.accumulate(a, src.to(dev), first=False, out=out)
    assert A.device_status() == A.FA_OK
    assert np.array_equal(a.cpu().numpy().view(np.uint32), want.view(np.uint32))
    assert torch.equal(out.cpu(), torch.from_numpy(want).to(torch.bfloat16))
    A.accumulate(a, src.to(dev), first=True)
    assert torch.equal(a.cpu(), src.float())
    out2 = torch.empty_like(out)
    A.accumulate(a, None, first=False, out=out2)                      # conversion only
    assert torch.equal(out2.cpu(), src) and torch.equal(a.cpu(), src.float())
    A.accumulate(a, None, first=True)                                 # zero
    assert not a.any()


def _problem(B, Hq, Hkv, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, h, N, D, generator=g).to(torch.bfloat16) for h in (Hq, Hkv, Hkv, Hq)]


def _virtual_ring(q, k, v, do, R, causal, scale):
    dev = _gpu()
    sh = lambda x: [cp.shard_sequence(x.to(dev), r, R) for r in range(R)]  # noqa: E731
    qs, ks, vs, dos = sh(q), sh(k), sh(v), sh(do)
    fw = cp.virtual_ring_fwd(qs, ks, vs, causal, scale)
    bw = cp.virtual_ring_bwd(qs, ks, vs, [f[0] for f in fw], dos, [f[1] for f in fw], causal, scale)
    assert A.device_status() == A.FA_OK, f"device status sites={A.timeout_sites():#x}"
    o = cp.unshard_sequence([f[0] for f in fw])
    lse = cp.unshard_sequence([f[1][..., None] for f in fw])[..., 0]
    grads = [cp.unshard_sequence([b[i] for b in bw]) for i in range(3)]
    return {n: _f64(t) for n, t in zip(("o", "lse", "dq", "dk", "dv"), [o, lse] + grads)}


CASES = [  # R, causal, B, Hq, Hkv, C, D
    (2, True, 1, 4, 2, 128, 128),
    (4, True, 1, 2, 2, 200, 64),      # chunks that are not a multiple of the 128-row tile
    (3, False, 2, 4, 1, 96, 128),
    (4, True, 1, 8, 8, 256, 128),
    (1, True, 1, 2, 1, 300, 128),     # one rank: the two chunks of the zigzag alone
]


@pytest.mark.parametrize("R,causal,B,Hq,Hkv,C,D", CASES)
def test_virtual_ring_matches_full_sequence(R, causal, B, Hq, Hkv, C, D):
    N = 2 * R * C
    q, k, v, do = _problem(B, Hq, Hkv, N, D, 1000 + R * 10 + D)
    scale = 1.0 / math.sqrt(D)
    g = _virtual_ring(q, k, v, do, R, causal, scale)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, scale, causal)
    dq_ref, dk_ref, dv_ref = oracle.attention_backward(q, k, v, do, scale, causal)
    assert np.abs(g["o"] - o_ref).max() <= O_TOL
    assert np.abs(g["lse"] - lse_ref).max() <= LSE_TOL
    for nm, ref in (("dq", dq_ref), ("dk", dk_ref), ("dv", dv_ref)):
        e = rel_fro(g[nm], ref)
        assert e <= G_TOL, f"{nm} rel Frobenius err {e}"


@pytest.mark.timeout(900)
def test_virtual_ring_long_sequence_sampled():
    """8 ranks' worth of a 16K-token GQA sequence (2048-row chunks), checked on
    sampled query and key rows of two K/V heads against the oracle."""
    R, B, Hq, Hkv, N, D = 4, 1, 8, 2, 16384, 128
    q, k, v, do = _problem(B, Hq, Hkv, N, D, 4242)
    scale = 1.0 / math.sqrt(D)
    g = _virtual_ring(q, k, v, do, R, True, scale)
    C = N // (2 * R)
    rows = np.array(sample_indices(N, 96, 9, must=(0, C - 1, C, 2 * C - 1, N // 2, N - C, N - 1)))
    for hkv in (0, 1):
        dq_s, dk_s, dv_s = oracle.attention_backward_sampled(q, k, v, do, scale, True, 0, hkv, rows, rows)
        G = Hq // Hkv
        for gi in range(G):
            h = hkv * G + gi
            o_r, lse_r = oracle.attention_forward_rows(q, k, v, scale, True, 0, h, rows)
            assert np.abs(g["o"][0, h, rows] - o_r).max() <= O_TOL
            assert np.abs(g["lse"][0, h, rows] - lse_r).max() <= LSE_TOL
            assert rel_fro(g["dq"][0, h, rows], dq_s[gi]) <= G_TOL
        assert rel_fro(g["dk"][0, hkv, rows], dk_s) <= G_TOL
        assert rel_fro(g["dv"][0, hkv, rows], dv_s) <= G_TOL
