"""float64 CPU arithmetic for the context-parallel schedule (tests only).

Plugs the oracle's per-pair forward, log-sum-exp merge and per-key-block
backward into tiled_attention_16_b200.context_parallel in place of the CUDA
kernels, so that the ring schedule, the zigzag layout and the exchange can be
checked on CPU (and over gloo) against the full-sequence oracle.
"""
import torch

import oracle


def _t(x):
    return torch.from_numpy(x)


class OracleOps:
    acc_dtype = torch.float64

    def empty_acc(self, shape, like):
        return torch.empty(shape, dtype=torch.float64, device=like.device)

    def fwd(self, q, k, v, causal_flag, scale):
        # a pair is either the causal diagonal (same positions) or entirely below it
        o, lse = oracle.attention_forward(q, k, v, scale, causal_flag)
        return _t(o), _t(lse)

    def bwd(self, q, k, v, o, do, lse, causal_flag, scale):
        dq, dk, dv = oracle.attention_backward_block(q, k, v, o, do, lse, scale, causal_flag, 0, 0)
        return _t(dq), _t(dk), _t(dv)

    def merge(self, o_acc, lse_acc, o_part, lse_part, first, out=None):
        if first:
            o_acc.copy_(o_part)
            lse_acc.copy_(lse_part)
        else:
            o, lse = oracle.merge_partials([o_acc, o_part], [lse_acc, lse_part])
            o_acc.copy_(_t(o))
            lse_acc.copy_(_t(lse))
        if out is not None:
            out.copy_(o_acc)

    def fwd_merge(self, q, k, v, causal_flag, scale, o_acc, lse_acc, first, out=None):
        o_p, lse_p = self.fwd(q, k, v, causal_flag, scale)
        self.merge(o_acc, lse_acc, o_p, lse_p, first, out)

    def bwd_prepare(self, o, do, lse, scale):
        # the oracle's block backward takes the full rows' output and LSE
        return (o, lse)

    def bwd_accumulate(self, q, k, v, do, prep, causal_flag, scale, dq_acc, dk_acc, dv_acc, first_dq, first_dkv):
        o, lse = prep
        dq, dk, dv = self.bwd(q, k, v, o, do, lse, causal_flag, scale)
        self.accumulate(dq_acc, dq, first_dq)
        self.accumulate(dk_acc, dk, first_dkv)
        self.accumulate(dv_acc, dv, first_dkv)

    def accumulate(self, acc, src, first, out=None):
        if first:
            acc.zero_()
        if src is not None:
            acc.add_(src)
        if out is not None:
            out.copy_(acc)
