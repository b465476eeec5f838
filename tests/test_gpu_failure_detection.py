"""Failure detection on the GPU, without a fault: a bounded wait that runs out.

fa_selftest_wait_timeout launches one CTA whose thread waits, with the same
bounded mbarrier wait every kernel of the library uses, on a barrier that
nothing completes.  After the wait limit (2 s) the wait must give up, record
its site in the device status word and raise the CTA abort flag; a second
waiter, started a quarter of the limit later, must leave through that flag
without recording its own site.  The host then reads FA_ERR_TIMEOUT with
exactly the first site, the word is cleared, and the context still computes
attention correctly.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    assert A.device_status(dev) == A.FA_OK          # nothing pending from earlier tests
    t0 = time.time()
    A.selftest_wait_timeout(site=5, site2=6)
    st = A.device_status(dev)                        # synchronises: the kernel ran about one wait limit
    waited = time.time() - t0
    assert st == A.FA_ERR_TIMEOUT
    assert A.timeout_sites() == 1 << 5               # the second waiter left through the abort flag
    assert 1.5 < waited < 60.0
    assert A.device_status(dev) == A.FA_OK           # the word was cleared
    # the context is still usable: a small forward against the oracle
    wl = Workload("after_timeout", B=1, Hq=2, Hkv=1, N=300, D=64, causal=True, seed=91)
    q, k, v, _ = make_inputs(wl)
    o, lse = A.fwd(q.to(dev), k.to(dev), v.to(dev), causal=True)
    assert A.device_status(dev) == A.FA_OK
    o_ref, lse_ref = oracle.attention_forward(q, k, v, wl.softmax_scale, True)
    assert np.abs(o.float().cpu().double().numpy() - o_ref).max() <= 2e-2
    assert np.abs(lse.double().cpu().numpy() - lse_ref).max() <= 1e-3
