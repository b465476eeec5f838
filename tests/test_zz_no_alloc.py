"""fa_bwd_noalloc: the backward entry point that allocates nothing.

Some callers cannot allocate device memory on the backward path: plugins whose
host runtime owns every device allocation, or latency-bound code where an
allocation is not acceptable.  fa_bwd_noalloc serves them with a fixed scratch
region the library reserves statically on each device.  This test calls it
through the C ABI twice in a row and checks each result against the regular
fa_bwd entry point (which takes a caller workspace) with the tolerance the
parity tests use.  The file is named to be collected last.
"""
import math

import numpy as np
import pytest
import torch

from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

G_TOL = 2e-2


def rel_fro(a, b):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * math.sqrt(b.size)))


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [(2, 8, 2, 1500, 128, True), (1, 4, 4, 333, 64, False)])
def test_noalloc_matches_workspace_backward_twice(B, Hq, Hkv, N, D, causal):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    wl = Workload("noalloc", B=B, Hq=Hq, Hkv=Hkv, N=N, D=D, causal=causal, seed=77)
    assert A.workspace_bytes(B, Hq, Hkv, N, D) <= A.NOALLOC_SCRATCH_BYTES
    q, k, v, do = (x.to(dev) for x in make_inputs(wl))
    o, lse = A.fwd(q, k, v, causal=causal)
    ref = A.bwd(q, k, v, o, do, lse, causal=causal)
    for call in range(2):
        got = A.bwd_noalloc(q, k, v, o, do, lse, causal=causal)
        assert A.device_status(dev) == A.FA_OK, f"call {call}: sites {A.timeout_sites():#x}"
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            e = rel_fro(g, r)
            assert e <= G_TOL, f"call {call}: {name} differs from fa_bwd, rel err {e}"


def test_noalloc_rejects_oversized_problem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    B, H, N, D = 1, 64, 81920, 64  # row statistics alone: 2 x 64 x 81920 x 4 B = 40 MiB
    assert A.workspace_bytes(B, H, H, N, D) > A.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(B, H, N, D, device=dev, dtype=torch.bfloat16)
    lse = torch.zeros(B, H, N, device=dev, dtype=torch.float32)
    with pytest.raises(A.FAError) as ei:
        A.bwd_noalloc(x, x, x, x, x, lse)
    assert ei.value.status == A.FA_ERR_TOO_LARGE
