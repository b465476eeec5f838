"""The kernels under CUDA-graph capture.

Launch-bound uses (small problems, one decode step per generated token) want
the launches captured once and replayed.  Every entry point enqueues only
kernels on the caller's stream and allocates nothing on the device, so a
forward + backward step and a decode call can be captured with
torch.cuda.graph and replayed.  In the deterministic backward mode each
replay must equal the eager result bit for bit, also after the inputs are
overwritten in place between replays; in the fused mode dQ is summed by fp32
reductions in varying order, so it is held to a tight relative error and
everything else to bitwise equality.
"""
import pytest
import torch

from tiled_attention_16_b200 import attention as A
from tiled_attention_16_b200.workloads import KvWorkload, Workload, make_inputs, make_kv_inputs

pytestmark = pytest.mark.gpu


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _rel(a, b):
    return float((a.float() - b.float()).norm() / b.float().norm().clamp_min(1e-6))


def _assert_replay(got_all, ref_all, fused):
    for i, (got, ref) in enumerate(zip(got_all, ref_all)):
        if fused and i == 2:   # dq
            assert _rel(got, ref) <= 2e-3
        else:
            assert torch.equal(got, ref)


@pytest.mark.parametrize("mode", ["deterministic", "fused"])
def test_forward_backward_step_replays(mode):
    dev = _gpu()
    with A.bwd_mode(mode):
        _step_replays(dev, mode == "fused")


def _step_replays(dev, fused):
    wl = Workload("graph", B=1, Hq=4, Hkv=2, N=1000, D=128, causal=True, seed=123)
    q, k, v, do = (x.to(dev) for x in make_inputs(wl))
    o, lse = torch.empty_like(q), torch.empty(1, 4, 1000, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(A.workspace_bytes(1, 4, 2, 1000, 128, True), device=dev, dtype=torch.uint8)

    def step():
        A.fwd(q, k, v, causal=True, out=o, lse=lse)
        A.bwd(q, k, v, o, do, lse, causal=True, dq=dq, dk=dk, dv=dv, workspace=ws)

    step()   # eager first: the library's one-time lookups happen outside capture
    torch.cuda.synchronize()
    eager = [t.clone() for t in (o, lse, dq, dk, dv)]
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream(dev).wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert A.device_status(dev) == A.FA_OK
    _assert_replay((o, lse, dq, dk, dv), eager, fused)
    # new inputs written in place: the replay computes on them
    q.copy_(torch.flip(q, dims=[2]))
    step()
    torch.cuda.synchronize()
    eager2 = [t.clone() for t in (o, lse, dq, dk, dv)]
    for t in (o, lse, dq, dk, dv):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert A.device_status(dev) == A.FA_OK
    _assert_replay((o, lse, dq, dk, dv), eager2, fused)
    assert not torch.equal(eager2[0], eager[0])


def test_decode_replays_bitwise():
    dev = _gpu()
    kw = KvWorkload("graph_kv", B=2, Hq=8, Hkv=2, Nq=1, Nk=5000, D=128, causal=True, seed=7)
    q, k, v = (x.to(dev) for x in make_kv_inputs(kw))
    o = torch.empty_like(q)
    lse = torch.empty(2, 8, 1, device=dev, dtype=torch.float32)
    ws = torch.empty(A.decode_workspace_bytes(2, 8, 2, 1, 5000, 128), device=dev, dtype=torch.uint8)

    def call():
        A.decode(q, k, v, causal=True, out=o, lse=lse, workspace=ws)

    call()
    torch.cuda.synchronize()
    ref_o, ref_l = o.clone(), lse.clone()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream(dev).wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    o.zero_()
    lse.zero_()
    for _ in range(5):
        g.replay()
    torch.cuda.synchronize()
    assert A.device_status(dev) == A.FA_OK
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)


def test_captured_forward_keeps_its_counter_slot():
    """A forward recorded into a CUDA graph takes a work-counter slot that no
    eager forward ever uses.  After more eager launches than the eager slot
    ring holds (so every eager slot has been reused), graph replays that run
    next to eager forwards on another stream still write every row, and both
    match their eager results bit for bit."""
    dev = _gpu()
    wl = Workload("graph_slot", B=2, Hq=8, Hkv=8, N=2048, D=128, causal=True, seed=31)
    q, k, v, _ = (x.to(dev) for x in make_inputs(wl))
    o_g = torch.empty_like(q)
    l_g = torch.empty(2, 8, 2048, device=dev, dtype=torch.float32)
    A.fwd(q, k, v, causal=True, out=o_g, lse=l_g)   # eager first: one-time lookups outside capture
    torch.cuda.synchronize()
    ref_o, ref_l = o_g.clone(), l_g.clone()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        A.fwd(q, k, v, causal=True, out=o_g, lse=l_g)
    torch.cuda.current_stream(dev).wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        A.fwd(q, k, v, causal=True, out=o_g, lse=l_g)
    torch.cuda.synchronize()
    # wrap the eager slot ring (1024 slots) with tiny forwards
    wt = Workload("tiny_slot", B=1, Hq=1, Hkv=1, N=128, D=64, causal=False, seed=32)
    tq, tk, tv, _ = (x.to(dev) for x in make_inputs(wt))
    for _ in range(1100):
        A.fwd(tq, tk, tv)
    torch.cuda.synchronize()
    # replays on one stream next to eager forwards of the same shape on another
    q2, k2, v2 = (torch.flip(x, dims=[2]).contiguous() for x in (q, k, v))
    ref2 = A.fwd(q2, k2, v2, causal=True)
    torch.cuda.synchronize()
    ref2 = tuple(t.clone() for t in ref2)
    side = torch.cuda.Stream(dev)
    outs = []
    for _ in range(6):
        o_g.zero_()
        l_g.zero_()
        torch.cuda.synchronize()
        g.replay()
        with torch.cuda.stream(side):
            for _ in range(4):
                outs.append(A.fwd(q2, k2, v2, causal=True))
        torch.cuda.synchronize()
        assert A.device_status(dev) == A.FA_OK
        assert torch.equal(o_g, ref_o) and torch.equal(l_g, ref_l)
    for o2, l2 in outs:
        assert torch.equal(o2, ref2[0]) and torch.equal(l2, ref2[1])
