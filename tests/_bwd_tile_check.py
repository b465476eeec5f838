"""Parity of the default (separate dQ pass) backward with the block of both
passes fixed by FA_BWD_TILE (m128: one CTA per 128 keys / query rows; m256: a
CTA pair per 256 keys / query rows with 256-row MMAs), run as a subprocess by test_gpu_parity.py because
the choice is read once per process.

Every case is compared with the fp64 oracle (relative Frobenius error of dQ,
dK, dV <= 2e-2); the list spans a pair whose second CTA has no keys, partial
key blocks in either CTA, the fully masked first query tile of the second
CTA, GQA/MQA groups and both masks.  Repeated calls must be bitwise equal.
Exits 0 when everything holds and the dK/dV and dQ kernels of the chosen block
ran, 1 otherwise.
"""
import math
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from tiled_attention_16_b200 import attention as A  # noqa: E402
from tiled_attention_16_b200.workloads import Workload, make_inputs  # noqa: E402

CASES = [  # B, Hq, Hkv, N, causal, sigma_qk
    (1, 2, 2, 1, True, 1.0), (1, 2, 1, 17, False, 1.0), (1, 2, 2, 128, True, 1.0), (1, 3, 3, 129, True, 1.0),
    (1, 4, 2, 200, True, 1.0), (2, 2, 2, 256, True, 1.0), (1, 4, 2, 257, False, 1.0), (1, 2, 2, 300, True, 3.0),
    (1, 8, 1, 384, True, 1.0), (1, 2, 2, 513, True, 1.0), (1, 4, 4, 640, False, 1.0), (1, 16, 2, 1000, True, 1.0),
    (2, 4, 2, 1500, True, 1.0),
]


def rel(g, r):
    g = g.float().cpu().double().numpy()
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-3 * math.sqrt(r.size)))


def main() -> int:
    tile = os.environ.get("FA_BWD_TILE", "")
    expect = {"m256": {"fa_bwd_dkdv_pair_kernel", "fa_bwd_dq_pair_kernel"},
              "m128": {"fa_bwd_dkdv_kernel", "fa_bwd_dq_kernel"}}[tile]
    dev = torch.device("cuda:0")
    A.set_bwd_mode("deterministic")   # the tile variants are those of the separate passes
    for (B, Hq, Hkv, N, causal, sqk) in CASES:
        wl = Workload("btile", B=B, Hq=Hq, Hkv=Hkv, N=N, D=128, causal=causal, seed=900 + N + Hq, sigma_qk=sqk)
        q, k, v, do = make_inputs(wl)
        sc = wl.softmax_scale
        qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
        o, lse = A.fwd(qd, kd, vd, causal=causal, scale=sc)
        A.profile_begin()
        g1 = A.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
        g2 = A.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
        ran = {name for name, (_, n) in A.profile_end().items() if n}
        if A.device_status(dev) != A.FA_OK or not expect <= ran:
            print(f"{tile}: bad status (sites {A.timeout_sites():#x}) or kernels {ran} for {wl}", flush=True)
            return 1
        if not all(torch.equal(a, b) for a, b in zip(g1, g2)):
            print(f"{tile}: repeated calls differ for {wl}", flush=True)
            return 1
        for name, g, r in zip(("dq", "dk", "dv"), g1, oracle.attention_backward(q, k, v, do, sc, causal)):
            e = rel(g, r)
            if e > 2e-2:
                print(f"{tile}: {name} rel err {e} for {wl}", flush=True)
                return 1
    print(f"{tile}: ok ({len(CASES)} shapes)", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
