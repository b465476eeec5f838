"""Parity of the backward in the dQ mode selected by FA_DQ_MODE (run as a
subprocess by test_gpu_parity.py; the mode is read once per process).

Exits 0 when every case matches the fp64 oracle within the parity tolerances
and the expected kernels ran, 1 otherwise.
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

CASES = [(1, 2, 2, 128, 64, False), (2, 3, 3, 17, 128, True), (1, 4, 2, 300, 128, True),
         (1, 8, 1, 384, 64, True), (1, 2, 2, 1, 128, True), (1, 16, 2, 256, 128, False)]


def main() -> int:
    mode = os.environ.get("FA_DQ_MODE", "auto")
    dev = torch.device("cuda:0")
    for (B, Hq, Hkv, N, D, causal) in CASES:
        wl = Workload("mode", B=B, Hq=Hq, Hkv=Hkv, N=N, D=D, causal=causal, seed=500 + N + D)
        q, k, v, do = make_inputs(wl)
        sc = wl.softmax_scale
        qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
        o, lse = A.fwd(qd, kd, vd, causal=causal, scale=sc)
        fused = mode in ("atomic", "fused") or (mode == "auto" and D == 128)   # auto: fused for D = 128
        expect = ({"fa_bwd_fused_kernel" if D == 128 else "fa_bwd_kernel", "fa_bwd_dq_convert"} if fused
                  else {"fa_bwd_dkdv_kernel", "fa_bwd_dq_kernel"})
        A.profile_begin()
        grads = A.bwd(qd, kd, vd, o, dod, lse, causal=causal, scale=sc)
        ran = {name for name, (_, n) in A.profile_end().items() if n}
        if A.device_status(dev) != A.FA_OK or not expect <= ran:
            print(f"{mode}: bad status or kernels {ran}", flush=True)
            return 1
        for name, g, r in zip(("dq", "dk", "dv"), grads, oracle.attention_backward(q, k, v, do, sc, causal)):
            g = g.float().cpu().double().numpy()
            e = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-3 * math.sqrt(r.size))
            if e > 2e-2:
                print(f"{mode}: {name} rel err {e} for {wl}", flush=True)
                return 1
    print(f"{mode}: ok", flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
