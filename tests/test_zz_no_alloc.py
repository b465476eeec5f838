"""fa_bwd_noalloc: the backward entry point that allocates nothing.

Some callers cannot allocate device memory on the backward path: plugins whose
host runtime owns every device allocation, or latency-bound code where an
allocation is not acceptable.  fa_bwd_noalloc serves them with a fixed scratch
region the library reserves statically on each device.  These tests call it
through the C ABI and check it:

  * twice in a row against the regular fa_bwd entry point (which takes a
    caller workspace) in its deterministic mode.  fa_bwd_noalloc always runs
    those passes, which have no floating-point reductions in global memory,
    so the two must agree bit for bit (unless FA_DQ_MODE forces the fused
    kernel on fa_bwd: then dQ, summed in varying order, is held to the parity
    tolerance instead);
  * once against the fp64 oracle at the parity tolerances;
  * after a call on a larger shape (ragged N, GQA, more rows of per-row
    statistics and a larger padded length) that leaves its contents in the
    shared scratch: the next, smaller call must still be exact.

The file is named to be collected last.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

G_TOL = 2e-2
FUSED = os.environ.get("FA_DQ_MODE") in ("atomic", "fused")   # the environment fixes fa_bwd's mode


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def rel_fro(a, b):
    a = a.float().cpu().double().numpy() if isinstance(a, torch.Tensor) else a
    b = b.float().cpu().double().numpy() if isinstance(b, torch.Tensor) else b
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-3 * math.sqrt(b.size)))


def assert_same(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        if FUSED and name == "dq":
            e = rel_fro(g, r)
            assert e <= G_TOL, f"{what}: {name} differs from fa_bwd, rel err {e}"
        else:
            assert torch.equal(g, r), f"{what}: {name} not bitwise equal to fa_bwd"


def inputs(dev, B, Hq, Hkv, N, D, causal, seed):
    wl = Workload("noalloc", B=B, Hq=Hq, Hkv=Hkv, N=N, D=D, causal=causal, seed=seed)
    with A.bwd_mode("deterministic"):   # the scratch fa_bwd_noalloc needs
        assert A.workspace_bytes(B, Hq, Hkv, N, D) <= A.NOALLOC_SCRATCH_BYTES
    cpu = make_inputs(wl)
    q, k, v, do = (x.to(dev) for x in cpu)
    o, lse = A.fwd(q, k, v, causal=causal)
    return cpu, (q, k, v, o, do, lse)


@pytest.mark.parametrize("B,Hq,Hkv,N,D,causal", [(2, 8, 2, 1500, 128, True), (1, 4, 4, 333, 64, False)])
def test_noalloc_matches_workspace_backward_twice(B, Hq, Hkv, N, D, causal):
    dev = _gpu()
    cpu, (q, k, v, o, do, lse) = inputs(dev, B, Hq, Hkv, N, D, causal, seed=77)
    with A.bwd_mode("deterministic"):
        ref = A.bwd(q, k, v, o, do, lse, causal=causal)
    for call in range(2):
        got = A.bwd_noalloc(q, k, v, o, do, lse, causal=causal)
        assert A.device_status(dev) == A.FA_OK, f"call {call}: sites {A.timeout_sites():#x}"
        assert_same(got, ref, f"call {call}")
    # and against the oracle (the exact gradients of the bf16 inputs)
    sc = 1.0 / math.sqrt(D)
    grads = oracle.attention_backward(cpu[0], cpu[1], cpu[2], cpu[3], sc, causal)
    for name, g, r in zip(("dq", "dk", "dv"), got, grads):
        e = rel_fro(g, r)
        assert e <= G_TOL, f"{name} vs oracle: rel err {e}"


def test_noalloc_after_larger_shape():
    """A larger call leaves its row statistics and counters in the shared
    scratch; a following smaller call (other padded length, other head count)
    must re-initialise what it reads and match fa_bwd exactly."""
    dev = _gpu()
    big = (2, 16, 4, 3001, 128, True)     # ragged N, GQA 4, Npad 3072
    small = (1, 3, 1, 257, 128, True)     # MQA, Npad 384, ragged last tile
    _, tb = inputs(dev, *big, seed=91)
    _, ts = inputs(dev, *small, seed=92)
    with A.bwd_mode("deterministic"):
        ref_small = A.bwd(*ts, causal=True)
        ref_big = A.bwd(*tb, causal=True)
    for rnd in range(2):
        got_big = A.bwd_noalloc(*tb, causal=True)
        got_small = A.bwd_noalloc(*ts, causal=True)
        assert A.device_status(dev) == A.FA_OK, f"round {rnd}: sites {A.timeout_sites():#x}"
        assert_same(got_big, ref_big, f"round {rnd}, larger shape")
        assert_same(got_small, ref_small, f"round {rnd}, smaller shape after the larger one")


def test_noalloc_rejects_oversized_problem():
    dev = _gpu()
    B, H, N, D = 1, 64, 81920, 64  # row statistics alone: 2 x 64 x 81920 x 4 B = 40 MiB
    with A.bwd_mode("deterministic"):
        assert A.workspace_bytes(B, H, H, N, D) > A.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(B, H, N, D, device=dev, dtype=torch.bfloat16)
    lse = torch.zeros(B, H, N, device=dev, dtype=torch.float32)
    with pytest.raises(A.FAError) as ei:
        A.bwd_noalloc(x, x, x, x, x, lse)
    assert ei.value.status == A.FA_ERR_TOO_LARGE
